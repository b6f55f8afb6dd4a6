#!/usr/bin/env python
"""Benchmark of the Fathom decode-step key scan on B200.

One step = the per-decode-step hot path over a resident bit-plane index:
plan (reverse water-filling) -> threshold pre-pass -> variable-depth
candidate scan -> radix top-k per query head -> union per KV head, for all
layer-head groups of the workload.  The index is built once (prefill,
``fathom_pack``) before timing; its build is timed separately and reported
under ``pack``.

Default workload: Qwen3-8B-shaped decode step at 1M tokens -- 36 layers x 8
KV heads = 288 groups, 128 channels, 4 query heads per group, 48 plane bits
per token, k = 512.  Keys, queries and sigma^2 are seeded synthetic data
(``long_context_decode_bit_b200.inputs``).  The 20.5 GB index is far larger
than L2, so no flush is needed between steps.

``--impl reference`` times the CPU oracle (test infrastructure) on the
host cores instead, on a bounded sample of the same workload.

Under torchrun every rank runs its own full workload (independent
sessions, weak scaling); only timing is reduced across ranks.
"""
from __future__ import annotations

import argparse
import dataclasses
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "keys scanned/s & scan GB/s vs HBM peak, 288 layer-heads @1M ctx, 48-bit"
FALLBACK_HBM_GBS = 6650.0


def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=("fathom", "reference"), default="fathom")
    ap.add_argument("--workload", default="qwen3-8b-step-288x1048576")
    ap.add_argument("--budget", type=int, default=48)
    ap.add_argument("--k", type=int, default=None)
    ap.add_argument("--no-sweep", action="store_true", help="skip the budget / per-layer sweep")
    ap.add_argument("--no-cpu", action="store_true", help="skip the CPU-oracle baseline")
    ap.add_argument("--cpu-groups", type=int, default=1, help="groups in the CPU-oracle sample")
    ap.add_argument("--host-resident", action="store_true",
                    help="index in page-locked host memory, read over the host link (multi-session case)")
    ap.add_argument("--sessions", type=int, default=3, help="sessions of the host-resident case")
    ap.add_argument("--case", choices=tuple(CASES), default=None,
                    help="one small timed case, for profiling a single kernel (see CASES)")
    ap.add_argument("--quiet", action="store_true")
    return ap.parse_args(argv)


# ----------------------------------------------------------------------------
# distributed plumbing (host logic; covered by tests with gloo on CPU)
# ----------------------------------------------------------------------------
def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", str(rank)))
    return rank, world, local


def rank_workload(w, rank: int):
    """Each rank scans its own independent sessions: same shapes, own seed."""
    return w if rank == 0 else dataclasses.replace(w, seed=w.seed + 7919 * rank)


def reduce_max(value: float, device=None) -> float:
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(device=None):
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        if device is not None and dist.get_backend() == "nccl":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


# ----------------------------------------------------------------------------
# clocks, peaks, profile-derived traffic
# ----------------------------------------------------------------------------
class ClockSampler:
    """nvidia-smi samples (every 50 ms) while the timed region runs."""
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.gpu_id = gpu_id
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.gpu_id, f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def _read(self):
        for ln in self.proc.stdout:
            self.lines.append(ln.strip())

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.thread.join(timeout=2)

    def summary(self):
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                smax = float(parts[1])
            except ValueError:
                continue
            for nm, v in zip(names, parts[4:8]):
                if v.lower().startswith("active"):
                    reasons.add(nm)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": smax, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": smax, "reasons": sorted(reasons),
                "samples": len(sm)}


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_HBM_GBS, "fallback"


def alu_roofline(fmas: int, ms: float, clocks: dict, props) -> dict:
    """The scan's binding roofline: its fp32 multiply-adds (G per key per
    active channel) against the FMA pipe, 128 lanes per SM per cycle at the
    SM clock sampled during the timed region."""
    mhz = clocks.get("sm_mhz") or clocks.get("sm_max_mhz") or 1965.0
    peak = props.multi_processor_count * 128 * mhz * 1e6 / 1e12
    achieved = fmas / (ms / 1e3) / 1e12
    return {"bound": "alu", "achieved": achieved, "peak": peak, "unit": "TFMA/s", "frac": achieved / peak,
            "what": "fp32 FMA pipe: SMs x 128 lanes x sampled SM clock; work = n x G x active channels",
            "fmas_per_launch": fmas}


def kernel_source_sha() -> str:
    h = hashlib.sha256()
    for name in ("scan.cu", "common.cuh", "ring.cuh"):
        with open(os.path.join(ROOT, "long_context_decode_bit_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def profiled_traffic(workload: str, budget: int):
    """DRAM bytes per launch of the filter scan from a committed ncu summary,
    if it was taken on the current kernel source; else None."""
    p = os.path.join(ROOT, "profiles", "scan_filter_traffic.json")
    try:
        with open(p) as f:
            d = json.load(f)
    except (OSError, ValueError):
        return None
    ent = d.get(f"{workload}@{budget}")
    if not ent or ent.get("kernel_sha") != kernel_source_sha():
        return None
    return float(ent["dram_bytes_per_launch"])


# ----------------------------------------------------------------------------
# GPU arm
# ----------------------------------------------------------------------------
def build_index(w, device, chunk: int = 8, log=print, rotated: bool = False):
    """Generate keys per chunk of groups and pack them at once (the raw keys
    of the full workload would not fit).  With ``rotated``, keys and
    queries are first expressed in each group's calibration eigenbasis.
    Returns planes, scales, sigma2, q and the pack timing of the second chunk."""
    import torch
    from long_context_decode_bit_b200 import basis, fathom, inputs
    nbs = fathom.nb_stride(w.n)
    planes = torch.zeros((w.H, w.D, 4, nbs), dtype=torch.int64, device=device)
    scales = torch.zeros((w.H, w.D, nbs), dtype=torch.int16, device=device)
    sigma2 = torch.empty((w.H, w.D), dtype=torch.float32, device=device)
    q = inputs.queries(w, 0, w.H, device=device).float().contiguous()
    pack_ms = None
    for h0 in range(0, w.H, chunk):
        h1 = min(w.H, h0 + chunk)
        keys = inputs.keys(w, h0, h1, device=device)
        U = None
        if rotated:
            # The basis and the rotated queries and calibration statistics are
            # small set-up work; the keys are rotated inside the pack kernel.
            U = basis.klt_basis(keys[:, :w.n_cal], q[h0:h1]).contiguous()
            q[h0:h1] = basis.rotate(q[h0:h1], U)
            sigma2[h0:h1] = inputs.calibration_sigma2(basis.rotate(keys[:, :w.n_cal], U), w.n_cal)
        else:
            sigma2[h0:h1] = inputs.calibration_sigma2(keys, w.n_cal)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        if rotated:
            fathom.pack_rotated(keys, U, planes=planes[h0:h1], scales=scales[h0:h1])
        else:
            fathom.pack(keys, planes=planes[h0:h1], scales=scales[h0:h1])
        e1.record()
        # Time the second chunk (the first launch of a kernel also loads it).
        if pack_ms is None and (h0 > 0 or h1 == w.H):
            torch.cuda.synchronize()
            pack_ms = (e0.elapsed_time(e1), h1 - h0, keys.numel() * keys.element_size())
        del keys
    torch.cuda.synchronize()
    ms, groups, kbytes = pack_ms
    out_bytes = groups * w.D * (4 * 8 + 2) * w.nb
    pack = {"ms_per_group": ms / groups, "keys_GBps": kbytes / ms / 1e6,
            "traffic_GBps": (kbytes + out_bytes) / ms / 1e6, "groups_timed": groups,
            "kernel": "pack_rotated_kernel (fused KLT rotation)" if rotated else "pack_kernel"}
    if rotated:   # D fused multiply-adds per coordinate per token
        pack["fma_T_per_s"] = groups * w.n * w.D * w.D / (ms / 1e3) / 1e12
    return planes, scales, sigma2, q, pack


def plan_bytes(step, w):
    """Algorithmic bytes of one filter scan: per group n*sum(t)/8 plane bytes,
    2 bytes per active channel per 64-token block, and the fp32 queries."""
    from long_context_decode_bit_b200 import accounting
    depth, _, n_active, _ = step.plan_out
    bits = depth.to("cpu").int().sum(dim=1).tolist()
    na = n_active.to("cpu").tolist()
    return accounting.step_scan_bytes(w.n, bits, na, w.G, w.D), bits, na


def time_steps(step_fn, steps, warmup, device, kernel_events=False):
    import torch
    for _ in range(warmup):
        step_fn(None)
    torch.cuda.synchronize(device)
    barrier(device)
    torch.cuda.synchronize(device)
    pairs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s0.record()
    for i in range(steps):
        step_fn(pairs[i])
    s1.record()
    torch.cuda.synchronize(device)
    total_ms = s0.elapsed_time(s1)
    kern_ms = [a.elapsed_time(b) for a, b in pairs] if kernel_events else []
    barrier(device)
    return total_ms, kern_ms


def run_gpu(args):
    import torch
    import torch.distributed as dist
    from long_context_decode_bit_b200 import fathom, inputs

    rank, world, local = dist_env()
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    log = (lambda *a: print(*a, file=sys.stderr, flush=True)) if (rank == 0 and not args.quiet) else (lambda *a: None)
    fathom.load()

    base = inputs.WORKLOADS[args.workload]
    if args.k is not None:
        base = dataclasses.replace(base, k=args.k)
    w = rank_workload(base, rank)
    B, k = args.budget, w.k
    t0 = time.time()
    planes, scales, sigma2, q, pack = build_index(w, device, log=log)
    log(f"[bench] index built in {time.time() - t0:.1f}s: {w.H} groups x {w.n} tokens, "
        f"{(planes.numel() * 8 + scales.numel() * 2) / 1e9:.2f} GB")

    step = fathom.Step(planes, scales, w.n, sigma2, w.G, k, budget=B)
    launches_per_step = 5   # plan, sample scan, tau, filter scan, top-k (the union runs inside it)

    def one(ev):
        step.run_plan(q)
        step.run_prepare(q)
        if ev is not None:
            ev[0].record()
        step.run_filter(q)
        if ev is not None:
            ev[1].record()
        step.run_topk()

    # Warm up once and make sure no group needs the dense rerun.
    one(None)
    torch.cuda.synchronize(device)
    fallback = step.repair(q)
    if fallback:
        log(f"[bench] {fallback} groups overflowed the candidate pass; their dense rerun is timed")

        def one(ev, _inner=one):  # noqa: F811
            _inner(ev)
            step.repair(q)

    alg_bytes, bits, na = plan_bytes(step, w)
    alg_fmas = w.n * w.G * sum(na)   # one fp32 multiply-add per (key, query head, active channel)
    props = torch.cuda.get_device_properties(device)
    gpu_id = f"GPU-{props.uuid}" if getattr(props, "uuid", None) else str(local)
    with ClockSampler(gpu_id) as clk:
        total_ms, filt_ms = time_steps(one, args.steps, args.warmup, device, kernel_events=True)
    clocks = clk.summary()
    idx, uni, cnt = step.topk_out
    bad_after = int((cnt < 0).sum().item())
    total_ms = reduce_max(total_ms, device)
    filt_mean = reduce_max(statistics.fmean(filt_ms), device)
    ms_per_step = total_ms / args.steps
    keys_per_step = world * w.H * w.n
    value = keys_per_step / (ms_per_step / 1e3)
    peak, peak_src = measured_peaks()
    achieved = alg_bytes / (filt_mean / 1e3) / 1e9
    traffic = profiled_traffic(base.name, B)

    # End to end through the public API: per step, queries H2D from pinned
    # host memory, the step, and its results D2H into pinned host memory.
    q_host = q.to("cpu").pin_memory()
    q_dev = torch.empty_like(q)
    res_host = [torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in step.topk_out]

    def e2e_step(_):
        q_dev.copy_(q_host, non_blocking=True)
        step.run_plan(q_dev)
        step.run_prepare(q_dev)
        step.run_filter(q_dev)
        step.run_topk()
        for hsrc, dev_t in zip(res_host, step.topk_out):
            hsrc.copy_(dev_t, non_blocking=True)
        torch.cuda.synchronize(device)
        if bool((res_host[2] < 0).any()):
            step.repair(q_dev)
            for hsrc, dev_t in zip(res_host, step.topk_out):
                hsrc.copy_(dev_t, non_blocking=True)
            torch.cuda.synchronize(device)

    e2e_ms, _ = time_steps(e2e_step, args.steps, max(3, args.warmup // 2), device)
    e2e_ms = reduce_max(e2e_ms, device) / args.steps
    h2d = q_host.numel() * q_host.element_size()
    d2h = sum(t.numel() * t.element_size() for t in res_host)

    sweep = None
    if not args.no_sweep and world == 1:   # the sweep is a single-GPU report; scaling runs time the step only
        sweep = run_sweep(w, planes, scales, sigma2, q, k, device, log)

    result = {
        "metric": METRIC, "value": value, "unit": "keys/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": {"workload": base.name, "layer_heads": w.H, "n": w.n, "head_dim": w.D, "gqa": w.G,
                   "budget_bits": B, "k": k, "key_dtype": "bf16", "basis": "raw",
                   "parallelism": "weak: independent sessions per GPU" if world > 1 else "single GPU",
                   "l2": "no flush: the 20 GB index is read once per step, far above the 126 MB L2"},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "traffic": traffic, "kernel": "scan_kernel<4> (FILTER)",
                     "peak_source": f"{peak_src} hbm_gbs (copy)"},
        "alu_roofline": alu_roofline(alg_fmas, filt_mean, clocks, props),
        "scan": {"ms": filt_mean, "GBps": achieved, "alg_bytes": alg_bytes,
                 "read_bits_per_token": alg_bytes * 8 / (w.H * w.n),
                 "plane_bits_mean": statistics.fmean(bits), "active_channels_mean": statistics.fmean(na),
                 "active_channels_range": [min(na), max(na)]},
        "e2e": {"value": keys_per_step / (e2e_ms / 1e3), "unit": "keys/s", "ms_per_step": e2e_ms,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": launches_per_step * args.steps + (3 * fallback * args.steps if fallback else 0),
        "clocks": clocks, "pack": pack, "fallback_groups": fallback, "overflow_after_timing": bad_after,
    }
    if sweep is not None:
        result["sweep"] = sweep
    if rank == 0 and not args.no_cpu:
        result["cpu_baseline"] = cpu_baseline(w, k, B, args.cpu_groups, device, log)
    if world > 1:
        dist.destroy_process_group()
    return result if rank == 0 else None


def h2d_bandwidth(device, nbytes=1 << 30, reps=10):
    """Best-of-10 pinned host -> device copy bandwidth (GB/s): the link roofline."""
    import torch
    src = torch.empty(nbytes, dtype=torch.uint8, pin_memory=True)
    dst = torch.empty(nbytes, dtype=torch.uint8, device=device)
    best = 0.0
    for _ in range(reps):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        dst.copy_(src, non_blocking=True)
        e1.record()
        torch.cuda.synchronize(device)
        best = max(best, nbytes / (e0.elapsed_time(e1) / 1e3) / 1e9)
    return best


def run_host_resident(args):
    """Multi-session decode step with every session's index in page-locked
    host memory, scanned zero-copy over the host link.  The pages' case is 16
    sessions of 256k..1M tokens (about 205 GB); the session count is scaled to
    the host's memory and reported."""
    import torch
    from long_context_decode_bit_b200 import fathom, inputs
    torch.cuda.set_device(0)
    device = torch.device("cuda", 0)
    log = (lambda *a: print(*a, file=sys.stderr, flush=True)) if not args.quiet else (lambda *a: None)
    fathom.load()
    lens = inputs.session_lengths(args.sessions, 262144, 1048576, seed=4242)
    sessions = []
    t0 = time.time()
    for si, n in enumerate(lens):
        w = inputs.Workload(f"session{si}", H=288, n=n, seed=500 + si)
        planes, scales, s2, q, _ = build_index(w, device, log=log)
        hp = torch.empty(planes.shape, dtype=planes.dtype, pin_memory=True)
        hs = torch.empty(scales.shape, dtype=scales.dtype, pin_memory=True)
        hp.copy_(planes)
        hs.copy_(scales)
        del planes, scales
        torch.cuda.empty_cache()
        sessions.append((w, hp, hs, s2, q))
    host_gb = sum(x[1].numel() * 8 + x[2].numel() * 2 for x in sessions) / 1e9
    log(f"[bench] {len(lens)} host-resident sessions {lens} ({host_gb:.1f} GB pinned) in {time.time() - t0:.0f}s")
    link = h2d_bandwidth(device)
    out = {}
    for name, kw in (("B48", dict(budget=48)), ("fixed136_r32", dict(fixed_r=32))):
        steps = [fathom.Step(hp, hs, w.n, s2, w.G, w.k, **kw) for (w, hp, hs, s2, q) in sessions]

        def one(ev):
            for st, (w, hp, hs, s2, q) in zip(steps, sessions):
                st.run(q, check_overflow=False)
        one(None)
        torch.cuda.synchronize(device)
        fb = sum(st.repair(q) for st, (w, _, _, _, q) in zip(steps, sessions))
        alg = sum(plan_bytes(st, w)[0] for st, (w, *_) in zip(steps, sessions))
        tot, _ = time_steps(one, args.steps, args.warmup, device)
        ms = tot / args.steps
        keys = sum(w.H * w.n for (w, *_) in sessions)
        out[name] = {"ms_per_step": ms, "keys_per_s": keys / (ms / 1e3), "alg_bytes": alg,
                     "link_GBps": alg / (ms / 1e3) / 1e9, "link_frac": alg / (ms / 1e3) / 1e9 / link,
                     "fallback_groups": fb}
        del steps
    return {"metric": "host-resident multi-session step: keys scanned/s and host-link GB/s vs measured H2D roofline",
            "value": out["B48"]["keys_per_s"], "unit": "keys/s", "n_gpus": 1, "steps": args.steps,
            "warmup": args.warmup, "higher_is_better": True, "dtype": "f32", "data": "synthetic",
            "config": {"workload": "host-resident sessions, Qwen3-8B shape (288 groups, D=128, G=4, k=512)",
                       "sessions": len(lens), "lengths": lens, "pinned_GB": host_gb,
                       "scaled_from": "16 sessions (about 205 GB) to fit the host's memory"},
            "link_roofline": {"h2d_GBps_best_of_10": link}, "budgets": out}


def run_sweep(w, planes, scales, sigma2, q, k, device, log):
    """Step time at other budgets, the fixed 136-bit scan on the same data,
    and the layer-sequential launch pattern (36 x 8 groups)."""
    import torch
    from long_context_decode_bit_b200 import fathom
    out = {}
    hbm_peak, _ = measured_peaks()
    fma_peak = torch.cuda.get_device_properties(device).multi_processor_count * 128 * 1965e6   # FMA lanes x max clock

    def fracs(moved_bytes, n, G, active, ms):
        """Filter scan's fraction of measured HBM bandwidth and of the fp32 FMA
        pipe (G multiply-adds per key per active channel, at the max SM clock)."""
        return {"hbm_frac": moved_bytes / (ms / 1e3) / 1e9 / hbm_peak,
                "fma_frac": n * G * sum(active) / (ms / 1e3) / fma_peak}
    variants = [(f"B{b}", dict(budget=b)) for b in (48, 68, 92, 136)] + [
        ("fixed136_r32", dict(fixed_r=32)),                        # 32 channels x 4 bits + scales
        ("sparq68_r16", dict(fixed_r=16)),                         # 16 channels x 4 bits + scales
        ("thumbnail_2bit", dict(fixed_r=w.D, fixed_bits=2))]       # 2 bits of every channel
    for name, kw in variants:
        st = fathom.Step(planes, scales, w.n, sigma2, w.G, k, **kw)

        def one(ev, st=st):
            st.run_plan(q)
            st.run_prepare(q)
            if ev is not None:
                ev[0].record()
            st.run_filter(q)
            if ev is not None:
                ev[1].record()
            st.run_topk()
        one(None)
        torch.cuda.synchronize(device)
        fb = st.repair(q)
        alg, bits, na = plan_bytes(st, w)
        tot, fk = time_steps(one, 5, 2, device, kernel_events=True)
        fm = statistics.fmean(fk)
        out[name] = {"ms_per_step": tot / 5, "scan_ms": fm, "scan_GBps": alg / (fm / 1e3) / 1e9,
                     "read_bits_per_token": alg * 8 / (w.H * w.n), "plane_bits_mean": statistics.fmean(bits),
                     "active_channels_mean": statistics.fmean(na), "fallback_groups": fb,
                     **fracs(alg, w.n, w.G, na, fm)}
        del st
    # The rotated-basis run on the Llama-3.1-8B shape (32 layers x 8 KV heads).
    from long_context_decode_bit_b200 import inputs as _inputs
    wl = _inputs.STEP_1M_LLAMA if w.n == _inputs.STEP_1M.n else dataclasses.replace(_inputs.STEP_1M_LLAMA, n=w.n)
    del_planes = None
    try:
        rp, rs, rs2, rq, rpack = build_index(wl, device, rotated=True)
        out["rotated_llama_pack"] = rpack
        for bname, bb in (("rotated_llama_B48", 48), ("rotated_llama_B136", 136)):
            st = fathom.Step(rp, rs, wl.n, rs2, wl.G, k, budget=bb)

            def one(ev, st=st):
                st.run_plan(rq)
                st.run_prepare(rq)
                if ev is not None:
                    ev[0].record()
                st.run_filter(rq)
                if ev is not None:
                    ev[1].record()
                st.run_topk()
            one(None)
            torch.cuda.synchronize(device)
            fb = st.repair(rq)
            alg, bits, na = plan_bytes(st, wl)
            tot, fk = time_steps(one, 5, 2, device, kernel_events=True)
            fm = statistics.fmean(fk)
            out[bname] = {"workload": wl.name, "ms_per_step": tot / 5, "scan_ms": fm,
                          "scan_GBps": alg / (fm / 1e3) / 1e9, "keys_per_s": wl.H * wl.n / (tot / 5 / 1e3),
                          "read_bits_per_token": alg * 8 / (wl.H * wl.n), "active_channels_mean": statistics.fmean(na),
                          "fallback_groups": fb, **fracs(alg, wl.n, wl.G, na, fm)}
            del st
        del rp, rs
        torch.cuda.empty_cache()
    except torch.cuda.OutOfMemoryError:
        out["rotated_llama"] = "skipped: not enough device memory"
    # Winner keys rebuilt from the planes for the union of the 48-bit step.
    st = fathom.Step(planes, scales, w.n, sigma2, w.G, k, budget=48)
    st.run(q)
    _, uni, cnt = st.topk_out
    rows_out = torch.empty((w.H, uni.shape[1], w.D), dtype=torch.float32, device=device)

    def rec(ev):
        fathom.dequant_rows(planes, scales, w.n, uni, cnt, out=rows_out)
    rec(None)
    tot, _ = time_steps(rec, 5, 2, device)
    nrows = int(cnt.clamp(min=0).sum().item())
    out["reconstruct_union_rows"] = {"ms": tot / 5, "rows": nrows, "rows_per_s": nrows / (tot / 5 / 1e3),
                                     "out_GBps": nrows * w.D * 4 / (tot / 5 / 1e3) / 1e9}
    # Per-layer budgets from the greedy split (mean 48 bits per group), on
    # the step's own queries and on an independent draw of calibration
    # queries, against the flat budget: step time and the relative expected
    # score error sum_l (sum_h sum_j w 4^-t / sum_h sum_j w) on the step's queries.
    from long_context_decode_bit_b200 import inputs as _inq
    nl = w.H // 8 if w.H % 8 == 0 else 1
    qf = q.float()
    wimp = sigma2 * (qf * qf).sum(1)

    def rel_err(budget):
        dp, _, _, _ = fathom.plan(sigma2, q, budget)
        e = (wimp.double() * torch.pow(4.0, -dp.double())).sum(1).view(nl, -1).sum(1)
        return float((e / wimp.double().sum(1).view(nl, -1).sum(1)).sum().item())
    q_cal = _inq.queries(dataclasses.replace(w, seed=w.seed + 1000), 0, w.H, device=device).float().contiguous()
    lb = {"layers": nl, "rel_error_flat": rel_err(48)}
    for tag, qc in (("in_sample", q), ("calibration_draw", q_cal)):
        bud = fathom.layer_budgets(sigma2, qc, nl, nl * 48)
        stl = fathom.Step(planes, scales, w.n, sigma2, w.G, k, budget=bud)

        def onel(ev, st=stl):
            st.run_plan(q)
            st.run_prepare(q)
            if ev is not None:
                ev[0].record()
            st.run_filter(q)
            if ev is not None:
                ev[1].record()
            st.run_topk()
        onel(None)
        torch.cuda.synchronize(device)
        fbl = stl.repair(q)
        tot, fk = time_steps(onel, 5, 2, device, kernel_events=True)
        bl = bud.view(nl, -1)[:, 0].tolist()
        lb[tag] = {"ms_per_step": tot / 5, "scan_ms": statistics.fmean(fk), "budget_min": min(bl),
                   "budget_max": max(bl), "rel_error": rel_err(bud), "fallback_groups": fbl}
        del stl
    out["per_layer_greedy_B48"] = lb
    # The fixed 136-bit scan over the nibble store (whole 4-bit codes): the
    # same bytes as the plane scan at depth 4, decoded from nibbles.
    nib = fathom.nibbles_from_planes(planes, w.n)
    stn = fathom.Step(planes, scales, w.n, sigma2, w.G, k, fixed_r=32, nibbles=nib)

    def onen(ev, st=stn):
        st.run_plan(q)
        st.run_prepare(q)
        if ev is not None:
            ev[0].record()
        st.run_filter(q)
        if ev is not None:
            ev[1].record()
        st.run_topk()
    onen(None)
    torch.cuda.synchronize(device)
    fbn = stn.repair(q)
    alg, bits, na = plan_bytes(stn, w)
    tot, fk = time_steps(onen, 5, 2, device, kernel_events=True)
    fm = statistics.fmean(fk)
    out["nibble136_r32"] = {"ms_per_step": tot / 5, "scan_ms": fm, "scan_GBps": alg / (fm / 1e3) / 1e9,
                            "read_bits_per_token": alg * 8 / (w.H * w.n), "fallback_groups": fbn,
                            **fracs(alg, w.n, w.G, na, fm)}
    del stn, nib
    torch.cuda.empty_cache()
    # The same scan over a token-major 4-bit copy (one D/2-byte row per token,
    # as a serving stack keeps a 4-bit K cache): whole rows move.
    from long_context_decode_bit_b200 import accounting as _acc
    tm = fathom.nibbles_tm_from_planes(planes, w.n)
    stt = fathom.Step(planes, scales, w.n, sigma2, w.G, k, fixed_r=32, nibbles=tm, token_major=True)

    def onet(ev, st=stt):
        st.run_plan(q)
        st.run_prepare(q)
        if ev is not None:
            ev[0].record()
        st.run_filter(q)
        if ev is not None:
            ev[1].record()
        st.run_topk()
    onet(None)
    torch.cuda.synchronize(device)
    fbt = stt.repair(q)
    na_t = stt.plan_out[2].to("cpu").tolist()
    alg_t = sum(_acc.token_major_scan_bytes(w.n, int(a), w.G, w.D) for a in na_t)
    useful = plan_bytes(stt, w)[0]
    tot, fk = time_steps(onet, 5, 2, device, kernel_events=True)
    fm = statistics.fmean(fk)
    out["nibble136_tm_r32"] = {"ms_per_step": tot / 5, "scan_ms": fm, "scan_GBps": alg_t / (fm / 1e3) / 1e9,
                               "moved_bits_per_token": alg_t * 8 / (w.H * w.n),
                               "useful_bits_per_token": useful * 8 / (w.H * w.n),
                               "store_bytes_per_token_per_kv_head": w.D // 2, "fallback_groups": fbt,
                               **fracs(alg_t, w.n, w.G, na_t, fm)}
    del stt, tm
    torch.cuda.empty_cache()
    # Attention of the step's query heads over their union rows, for the
    # first layer's 8 groups (their full-precision K/V cache regenerated).
    from long_context_decode_bit_b200 import inputs as _inp
    la = min(8, w.H)
    kc = _inp.keys(w, 0, la, device=device)
    vc = _inp.values(w, 0, la, device=device)
    uni8, cnt8 = uni[:la].contiguous(), cnt[:la].contiguous()
    q8 = q[:la].float().contiguous()
    att_out = torch.empty((la, w.G, w.D), dtype=torch.float32, device=device)
    att_ws = torch.empty(fathom.union_attention_workspace_bytes(la, w.G, w.D, uni8.shape[1]), dtype=torch.uint8,
                         device=device)

    def att(ev):
        fathom.union_attention(kc, vc, q8, uni8, cnt8, out=att_out, workspace=att_ws)
    att(None)
    tot, _ = time_steps(att, 5, 2, device)
    arows = int(cnt8.clamp(min=0).sum().item())
    out["union_attention_one_layer"] = {"groups": la, "ms": tot / 5, "rows": arows,
                                        "kv_bytes": arows * 2 * w.D * kc.element_size(),
                                        "kv_GBps": arows * 2 * w.D * kc.element_size() / (tot / 5 / 1e3) / 1e9}
    # The same kernel across a whole step's 288 groups: a 131,072-key K/V
    # cache per group and 2,048 scattered union rows each (random, sorted).
    aw = dataclasses.replace(w, name="attention-288x131072", n=131072, seed=w.seed + 7)
    try:
        kc2 = _inp.keys(aw, 0, aw.H, device=device)
        vc2 = _inp.values(aw, 0, aw.H, device=device)
        gen = torch.Generator(device=device)
        gen.manual_seed(97)
        M2 = w.G * k
        uni2 = torch.sort(torch.randperm(aw.n, generator=gen, device=device)[:M2].repeat(aw.H, 1), dim=1)[0]
        uni2 = uni2.to(torch.int32).contiguous()
        cnt2 = torch.full((aw.H,), M2, dtype=torch.int32, device=device)
        out2 = torch.empty((aw.H, w.G, w.D), dtype=torch.float32, device=device)
        ws2 = torch.empty(fathom.union_attention_workspace_bytes(aw.H, w.G, w.D, M2), dtype=torch.uint8, device=device)

        q2 = q.float().contiguous()

        def att2(ev):
            fathom.union_attention(kc2, vc2, q2, uni2, cnt2, out=out2, workspace=ws2)
        att2(None)
        tot, _ = time_steps(att2, 5, 2, device)
        nb2 = aw.H * M2 * 2 * w.D * kc2.element_size()
        out["union_attention_288_groups"] = {"groups": aw.H, "n": aw.n, "rows_per_group": M2, "ms": tot / 5,
                                             "kv_bytes": nb2, "kv_GBps": nb2 / (tot / 5 / 1e3) / 1e9}
        del kc2, vc2, uni2, cnt2, out2, ws2, q2
    except torch.cuda.OutOfMemoryError:
        out["union_attention_288_groups"] = "skipped: not enough device memory"
    del st, rows_out, kc, vc, att_out, att_ws
    # Session calibration from the session's own keys: one layer's 8 KV heads
    # and one KV head at n = 100,000, with and without the covariance.
    from long_context_decode_bit_b200 import inputs as _inputs
    cw = dataclasses.replace(_inputs.STEP_1M, name="calibration-8x100000", H=8, n=100_000, seed=21)
    ck = _inputs.keys(cw, 0, cw.H, device=device)
    cws = torch.empty(fathom.calibrate_workspace_bytes(cw.H, cw.D, True), dtype=torch.uint8, device=device)
    cal = {}
    for label, kk, cov in (("layer_8_heads_cov", ck, True), ("layer_8_heads_sigma2", ck, False),
                           ("one_head_cov", ck[:1], True)):
        def calf(ev, kk=kk, cov=cov):
            fathom.calibrate(kk, with_cov=cov, workspace=cws)
        calf(None)
        tot, _ = time_steps(calf, 5, 2, device)
        cal[label] = {"ms": tot / 5, "heads": kk.shape[0], "n": cw.n}
    out["calibrate_100k"] = cal
    del ck, cws
    layers = w.H // 8 if w.H % 8 == 0 else 1
    per = w.H // layers
    steps = [fathom.Step(planes[l * per:(l + 1) * per], scales[l * per:(l + 1) * per], w.n,
                         sigma2[l * per:(l + 1) * per], w.G, k, budget=48) for l in range(layers)]
    qs = [q[l * per:(l + 1) * per] for l in range(layers)]

    def seq(ev):
        for st, ql in zip(steps, qs):
            st.run(ql, check_overflow=False)
    seq(None)
    tot, _ = time_steps(seq, 5, 2, device)
    # The same launches replayed from a CUDA graph (no host issue cost).
    side = torch.cuda.Stream(device)
    side.wait_stream(torch.cuda.current_stream(device))
    with torch.cuda.stream(side):
        seq(None)
    torch.cuda.current_stream(device).wait_stream(side)
    torch.cuda.synchronize(device)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        seq(None)
    tg, _ = time_steps(lambda ev: graph.replay(), 5, 2, device)
    del graph
    out["per_layer_B48"] = {"layers": layers, "groups_per_layer": per, "ms_per_step": tot / 5,
                            "ms_per_step_graph": tg / 5, "launches_per_layer": 5}
    del steps
    out["host_resident_1M"] = host_resident_entry(w, planes, scales, sigma2, q, k, device, log)
    return out


def host_resident_entry(w, planes, scales, sigma2, q, k, device, log):
    """One session of the step's index (288 groups x 2^20 tokens, about 20 GB)
    in page-locked host memory, scanned zero-copy over the host link at B = 48
    and B = 136; bytes read per step against the measured H2D bandwidth
    (best of 10), with the clocks of the timed region."""
    import torch
    from long_context_decode_bit_b200 import fathom
    t0 = time.time()
    hp = torch.empty(planes.shape, dtype=planes.dtype, pin_memory=True)
    hs = torch.empty(scales.shape, dtype=scales.dtype, pin_memory=True)
    hp.copy_(planes)
    hs.copy_(scales)
    pinned_gb = (hp.numel() * 8 + hs.numel() * 2) / 1e9
    log(f"[bench] host-resident session: {pinned_gb:.1f} GB pinned in {time.time() - t0:.0f}s")
    link = h2d_bandwidth(device)
    props = torch.cuda.get_device_properties(device)
    gpu_id = f"GPU-{props.uuid}" if getattr(props, "uuid", None) else str(device.index or 0)
    out = {"workload": w.name, "pinned_GB": pinned_gb, "h2d_GBps_best_of_10": link}
    for bname, bb in (("B48", 48), ("B136", 136)):
        st = fathom.Step(hp, hs, w.n, sigma2, w.G, k, budget=bb)

        def one(ev, st=st):
            st.run(q, check_overflow=False)
        one(None)
        torch.cuda.synchronize(device)
        fb = st.repair(q)
        alg = plan_bytes(st, w)[0]
        with ClockSampler(gpu_id) as clk:
            tot, _ = time_steps(one, 6, 1, device)
        ms = tot / 6
        out[bname] = {"ms_per_step": ms, "keys_per_s": w.H * w.n / (ms / 1e3), "alg_bytes": alg,
                      "read_bits_per_token": alg * 8 / (w.H * w.n), "link_GBps": alg / (ms / 1e3) / 1e9,
                      "link_frac": alg / (ms / 1e3) / 1e9 / link, "fallback_groups": fb, "clocks": clk.summary()}
        del st
    del hp, hs
    return out


# ----------------------------------------------------------------------------
# CPU oracle (baseline leg and reference arm)
# ----------------------------------------------------------------------------
def _oracle_sample(w, groups: int, device):
    import numpy as np
    import torch
    import oracle
    from long_context_decode_bit_b200 import inputs
    k = inputs.keys(w, 0, groups, device=device)
    s2 = inputs.calibration_sigma2(k, w.n_cal).cpu().numpy()
    qn = inputs.queries(w, 0, groups, device=device).float().cpu().numpy()
    kn = k.contiguous().view(torch.int16).cpu().numpy().view(np.uint16) if k.dtype == torch.bfloat16 \
        else k.cpu().numpy()
    del k
    planes, scales = oracle.pack(kn)
    return planes, scales, s2, qn


def _oracle_step(planes, scales, s2, qn, n, B, k):
    import oracle
    depth = oracle.plan(s2, qn, B)[0]
    sc = oracle.scan(planes, scales, depth, qn, n, with_l1=False)
    oracle.topk(sc, k)


def _cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for ln in f:
                if ln.startswith("model name"):
                    return ln.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def _oracle_group_worker(args):
    """One process: oracle pack (untimed), then plan + scan + top-k of one group (timed)."""
    wname, seed, h, B, k = args
    import numpy as np
    import torch
    import oracle
    from long_context_decode_bit_b200 import inputs
    torch.set_num_threads(1)
    w = dataclasses.replace(inputs.WORKLOADS[wname], seed=seed)
    kk = inputs.keys(w, h, h + 1)
    s2 = inputs.calibration_sigma2(kk, w.n_cal).numpy()
    qn = inputs.queries(w, h, h + 1).float().numpy()
    kn = kk.contiguous().view(torch.int16).numpy().view(np.uint16) if kk.dtype == torch.bfloat16 else kk.numpy()
    planes, scales = oracle.pack(kn)
    t = time.perf_counter()
    _oracle_step(planes, scales, s2, qn, w.n, B, k)
    return time.perf_counter() - t


def cpu_baseline(w, k, B, groups, device, log):
    """The oracle on the host cores: one group on one core, then one group
    per core on every core at once (independent groups, separate processes)."""
    import multiprocessing as mpr
    planes, scales, s2, qn = _oracle_sample(w, groups, device)
    t = time.perf_counter()
    _oracle_step(planes, scales, s2, qn, w.n, B, k)
    dt = time.perf_counter() - t
    one_core = groups * w.n / dt
    cores = os.cpu_count() or 1
    all_cores = None
    try:
        ctx = mpr.get_context("spawn")
        jobs = [(w.name, w.seed, h, B, k) for h in range(min(cores, w.H))]
        t = time.perf_counter()
        with ctx.Pool(len(jobs)) as pool:
            times = pool.map(_oracle_group_worker, jobs)
        wall = time.perf_counter() - t
        all_cores = len(jobs) * w.n / max(times)   # slowest process bounds the parallel rate
        log(f"[bench] CPU oracle: 1 core {one_core / 1e6:.2f} M keys/s; {len(jobs)} cores "
            f"{all_cores / 1e6:.2f} M keys/s (wall incl. set-up {wall:.0f}s)")
    except Exception as e:   # a pool failure must not cost the GPU measurement
        log(f"[bench] all-core oracle run failed: {e}")
    use_all = all_cores is not None
    return {"value": all_cores if use_all else one_core, "unit": "keys/s",
            "cores": min(cores, w.H) if use_all else 1, "kind": "oracle",
            "single_core_value": one_core, "cpu_model": _cpu_model(), "nproc": cores,
            "sample": (f"plan + fp64 scan + full-sort top-k + union of whole groups at full length n={w.n} "
                       f"(keys packed by the oracle outside the timed region): one group per process on "
                       f"{min(cores, w.H)} processes at once, rate bounded by the slowest; single-core: "
                       f"{groups} group(s) on one core")}


def reference_keys(n: int, steps: int, warmup: int, groups: int, budget_s: float = 120.0,
                   keys_per_s: float = 0.6e6) -> int:
    """Keys per group of one reference-arm step: all n, or a prefix (whole
    2,048-key tiles, at least 8 of them) small enough that steps + warmup
    steps of the single-core oracle (about 0.6 M keys/s) take about budget_s."""
    n_s = int(budget_s * keys_per_s / max(1, steps + warmup) / max(1, groups)) // 2048 * 2048
    return max(min(n, n_s), min(n, 8 * 2048))


def run_reference(args):
    import torch
    rank, world, _ = dist_env()
    if rank != 0:
        return None
    from long_context_decode_bit_b200 import inputs
    base = inputs.WORKLOADS[args.workload]
    if args.k is not None:
        base = dataclasses.replace(base, k=args.k)
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    groups = max(1, args.cpu_groups)
    n_s = reference_keys(base.n, args.steps, args.warmup, groups)
    wl = dataclasses.replace(base, n=n_s) if n_s < base.n else base
    planes, scales, s2, qn = _oracle_sample(wl, groups, dev)
    for _ in range(args.warmup):
        _oracle_step(planes, scales, s2, qn, wl.n, args.budget, base.k)
    t = time.perf_counter()
    for _ in range(args.steps):
        _oracle_step(planes, scales, s2, qn, wl.n, args.budget, base.k)
    dt = (time.perf_counter() - t) / args.steps
    value = groups * wl.n / dt
    sample = (f"each step: {groups} of {base.H} groups, their first {wl.n} of n={base.n} keys (plan + fp64 scan + "
              f"full-sort top-k + union), single-threaded C oracle")
    return {"impl": "reference", "metric": METRIC, "value": value, "unit": "keys/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": base.name, "layer_heads": base.H, "n": base.n, "head_dim": base.D,
                       "gqa": base.G, "budget_bits": args.budget, "k": base.k},
            "cpu_baseline": {"value": value, "unit": "keys/s", "cores": 1, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "keys/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


# ----------------------------------------------------------------------------
# Small single-kernel cases (profiling targets; a few GB on the device)
# ----------------------------------------------------------------------------
def _case_layer(args, dev):
    """One layer of the step: 8 groups x 2^20 keys, B = 48 (the chain the
    layer-sequential step launches 36 times)."""
    from long_context_decode_bit_b200 import fathom, inputs
    w = dataclasses.replace(inputs.STEP_1M, H=8)
    planes, scales, s2, q, _ = build_index(w, dev, log=lambda *a: None)
    st = fathom.Step(planes, scales, w.n, s2, w.G, w.k, budget=48)
    return w, (lambda ev: st.run(q, check_overflow=False))


def _case_rows(args, dev):
    """The union's winner rows rebuilt from the planes, 288 groups x 131,072 keys."""
    import torch
    from long_context_decode_bit_b200 import fathom, inputs
    w = inputs.STEP_128K
    planes, scales, s2, q, _ = build_index(w, dev, log=lambda *a: None)
    st = fathom.Step(planes, scales, w.n, s2, w.G, w.k, budget=48)
    st.run(q)
    _, uni, cnt = st.topk_out
    out = torch.empty((w.H, uni.shape[1], w.D), dtype=torch.float32, device=dev)
    return w, (lambda ev: fathom.dequant_rows(planes, scales, w.n, uni, cnt, out=out))


def _case_attention(args, dev):
    """Attention over 2,048 scattered union rows per group, 32 groups of a
    131,072-key bf16 K/V cache."""
    import torch
    from long_context_decode_bit_b200 import fathom, inputs
    w = dataclasses.replace(inputs.STEP_1M, name="attention-32x131072", H=32, n=131072, seed=inputs.STEP_1M.seed + 7)
    kc, vc = inputs.keys(w, 0, w.H, device=dev), inputs.values(w, 0, w.H, device=dev)
    q = inputs.queries(w, 0, w.H, device=dev).float().contiguous()
    gen = torch.Generator(device=dev)
    gen.manual_seed(97)
    M = w.G * w.k
    uni = torch.sort(torch.randperm(w.n, generator=gen, device=dev)[:M].repeat(w.H, 1), dim=1)[0].to(torch.int32)
    cnt = torch.full((w.H,), M, dtype=torch.int32, device=dev)
    out = torch.empty((w.H, w.G, w.D), dtype=torch.float32, device=dev)
    ws = torch.empty(fathom.union_attention_workspace_bytes(w.H, w.G, w.D, M), dtype=torch.uint8, device=dev)
    return w, (lambda ev: fathom.union_attention(kc, vc, q, uni.contiguous(), cnt, out=out, workspace=ws))


def _case_token_major(args, dev):
    """The fixed 136-bit step over the token-major 4-bit copy, 16 groups x 2^20 keys."""
    from long_context_decode_bit_b200 import fathom, inputs
    w = dataclasses.replace(inputs.STEP_1M, H=16)
    planes, scales, s2, q, _ = build_index(w, dev, log=lambda *a: None)
    tm = fathom.nibbles_tm_from_planes(planes, w.n)
    st = fathom.Step(planes, scales, w.n, s2, w.G, w.k, fixed_r=32, nibbles=tm, token_major=True)
    return w, (lambda ev: st.run(q, check_overflow=False))


def _case_pack_rotated(args, dev):
    """Keys rotated inside the pack kernel: 8 Llama-shaped groups x 2^20 bf16 keys."""
    import torch
    from long_context_decode_bit_b200 import basis, fathom, inputs
    w = dataclasses.replace(inputs.STEP_1M_LLAMA, H=8)
    keys = inputs.keys(w, 0, w.H, device=dev)
    q = inputs.queries(w, 0, w.H, device=dev).float().contiguous()
    U = basis.klt_basis(keys[:, :w.n_cal], q).contiguous()
    nbs = fathom.nb_stride(w.n)
    planes = torch.zeros((w.H, w.D, 4, nbs), dtype=torch.int64, device=dev)
    scales = torch.zeros((w.H, w.D, nbs), dtype=torch.int16, device=dev)
    return w, (lambda ev: fathom.pack_rotated(keys, U, planes=planes, scales=scales))


CASES = {"pack-rotated-8x1048576": _case_pack_rotated, "layer-8x1048576": _case_layer, "rows-288x131072": _case_rows, "attention-32x131072": _case_attention,
         "token-major-16x1048576": _case_token_major}


def run_case(args):
    import torch
    from long_context_decode_bit_b200 import fathom
    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    fathom.load()
    w, fn = CASES[args.case](args, dev)
    fn(None)
    torch.cuda.synchronize(dev)
    tot, _ = time_steps(fn, args.steps, args.warmup, dev)
    return {"case": args.case, "workload": w.name, "steps": args.steps, "warmup": args.warmup,
            "ms_per_call": tot / args.steps}


def main(argv=None):
    args = parse_args(argv)
    if args.case is not None:
        res = run_case(args)
    elif args.impl == "reference":
        res = run_reference(args)
    elif args.host_resident:
        res = run_host_resident(args)
    else:
        res = run_gpu(args)
    if res is not None:
        print(json.dumps(res), flush=True)


if __name__ == "__main__":
    main()
